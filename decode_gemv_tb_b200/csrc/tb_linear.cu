// tb_linear.cu -- y = W x (and Y = X W^T for M <= 16) straight from the
// packed 2- and 3-bit codewords.
//
// ThinkBit page "ThinkBit은 2비트 양자화에서 추론 능력 보존을 추론 평가로
// 검증한다" (onedev.kr/papers/1416): section 무엇인가 -- every decoded token
// reads every weight, so decode is bound by memory bandwidth; section
// 어떻게 동작하나 -- w = c * s, one bf16 scale per 128 weights, dequant is one
// multiply; section 전제와 한계 -- no kernel read the 2/3-bit codes directly,
// which is why checkpoints ship in 4-bit containers.
//
// The arithmetic per output row n and 128-group g is
//     y[n] += s[n][g] * (sum_k u[n][k] x[k]  -  offset * sum_k x[k])
// with u = c + offset the stored code (offset 2 or 4), so the codes never
// need to be turned into signed values; the second sum does not depend on
// the row and is computed once per call.
//
// Decode without arithmetic.  A bf16 bit pattern P < 256 (exponent field 0
// or 1) has the value P * 2^-133 exactly.  Masking one 2-bit field at bit
// position p of each 16-bit half of a packed word therefore yields a bf16x2
// register holding u * 2^(p-133) for two codes: one LOP3 per code pair, no
// conversion, no magic-number subtraction.  The factor 2^(133-p) is folded
// into the activations: a small preparation kernel writes
//     xs[k] = x[k] * 2^(133 - S_g - p(k))          (exact: powers of two)
// where S_g = exponent(max |x| of group g) + 7 keeps xs inside the bf16
// range, plus per group (offset * sum x, 2^S_g).  The tensor pipe then
// computes sum u * x * 2^-S_g exactly product by product, accumulating in
// fp32 (mma.sync m16n8k16 bf16, the multiply-accumulate off the ALU and FMA
// pipes, which the decode needs: at 2.125 bits/weight the SM has about 0.7
// integer-pipe operations per weight at full HBM speed).
//
// Work split: a CTA of 8 warps owns 8/S tiles of 16 rows; the S warps of a
// tile split K by contiguous 128-groups and reduce through shared memory in
// a fixed order (deterministic, no atomics, no scratch beyond the prepared
// activations).  Each warp streams its rows' packed codes into a private
// shared-memory ring with L1-bypassing cp.async copies, kStages - 1 groups
// ahead, so no registers are held by loads in flight.  The main kernel is a
// programmatic dependent of the preparation kernel: it starts its weight
// copies before waiting for the prepared activations.
#include "tb_device.cuh"
#include "tb_internal.h"
#include "tb_partition.h"

#include <algorithm>

namespace tb {
namespace {

constexpr int kWarps = 8;
constexpr int kThreads = kWarps * 32;

// ---- decode tables ---------------------------------------------------------
// A decoded register holds the stored codes u of two codes as
// bf16 u * 2^(p - 133): p is the field's bit position inside its 16-bit half
// after masking.  The preparation kernel multiplies each activation by
// 2^(133 - S - p) of the field its code lands in, and stores the activations
// in the order the MMAs consume them.
//
// 2-bit word (16 codes k = 0..15, field m = codes 2m, 2m+1 at bits 2m and
// 16+2m): fields 0..3 masked in place (p = 2m), fields 4..7 after >> 8
// (p = 2m - 8).  MMA r of a word takes fields 2r, 2r+1 = codes 4r .. 4r+3,
// natural order.
__device__ __forceinline__ int pos_int2(int m) { return 2 * (m & 3); }

// 3-bit block (32 codes, field m = codes 2m, 2m+1 = bit m / 16+m of each
// plane).  Field positions after the decode below, and the two fields each
// of the eight MMAs takes (A-operand k-slots 0-1 and 8-9 hold the first
// field, 2-3 and 10-11... i.e. register a0/a1 = first field, a2/a3 = second).
__constant__ int8_t kPosInt3[16] = {0, 1, 2, 3, 4, 5, 0, 1, 2, 3, 4, 5, 0, 1, 0, 1};
__constant__ int8_t kMmaFieldInt3[8][2] = {{0, 1}, {3, 4}, {6, 7}, {9, 10}, {12, 13}, {2, 5}, {8, 11}, {14, 15}};

__device__ __forceinline__ uint32_t shr_fma(uint32_t x, int k) { return __umulhi(x, 1u << (32 - k)); }

// masks with a bit at first + 3i + shift (i < count) in both halves
constexpr uint32_t bits_at(int first, int count, int shift) {
    uint32_t m = 0;
    for (int i = 0; i < count; ++i) m |= (1u << (first + 3 * i + shift)) | (1u << (16 + first + 3 * i + shift));
    return m;
}

// d = A B (first MMA of a group: C is the constant zero, no re-zeroing of d)
__device__ __forceinline__ void mma16816_z(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                           uint32_t b0, uint32_t b1) {
    asm volatile(
        "{\n .reg .f32 z;\n mov.f32 z, 0f00000000;\n"
        " mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {z,z,z,z};\n}"
        : "=f"(d[0]), "=f"(d[1]), "=f"(d[2]), "=f"(d[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

__device__ __forceinline__ void mma16816(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                         uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%0,%1,%2,%3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// ---- cp.async (global -> shared, L1 bypass) ---------------------------------------
__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(dst), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_wait() {
    asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}
__device__ __forceinline__ uint32_t smem_u32(const void* p) { return (uint32_t)__cvta_generic_to_shared(p); }

// ---------------------------------------------------------------------------
// Preparation: one warp per (item, activation row m, group g).
__global__ void __launch_bounds__(kThreads) k_prep(const __grid_constant__ Launch L, int total_warps) {
    pdl_trigger();  // the main kernel may start streaming weights now
    const int wi = blockIdx.x * kWarps + (threadIdx.x >> 5), lane = threadIdx.x & 31;
    if (L.zero) {  // stream-K tile counters (the previous call may still use them: after the wait)
        pdl_wait();
        for (int i = blockIdx.x * kThreads + threadIdx.x; i < L.n_zero; i += gridDim.x * kThreads) L.zero[i] = 0;
    }
    if (wi >= total_warps) return;
    int ii = 0;
    for (int i = 1; i < L.n_items; ++i)
        if (wi >= L.it[i].prep_begin) ii = i;
    const Item& I = L.it[ii];
    const int64_t K = I.K;
    const int M = I.M, grid = I.grid;
    const int64_t wl = wi - I.prep_begin;
    const int64_t grp = wl / M;
    const int m = (int)(wl - grp * M);
    pdl_wait();  // x may be written by the previous kernel in the stream
    const uint16_t* xg = I.X + m * I.ldx + grp * kGroup;
    // group statistics over the natural order: lane holds x[4 lane .. 4 lane + 3]
    const uint2 raw = __ldg(reinterpret_cast<const uint2*>(xg + 4 * lane));
    const uint32_t hv[4] = {raw.x & 0xFFFFu, raw.x >> 16, raw.y & 0xFFFFu, raw.y >> 16};
    int e = 0;
    float sum = 0.f;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        e = max(e, (int)((hv[j] >> 7) & 0xFFu));
        sum += bf16_bits_to_float(hv[j]);
    }
#pragma unroll
    for (int o = 16; o; o >>= 1) {
        e = max(e, __shfl_xor_sync(0xffffffffu, e, o));
        sum += __shfl_xor_sync(0xffffffffu, sum, o);
    }
    // S = exponent of max|x| + 7 (a zero / subnormal group counts as 2^-126)
    const int S = min(max(e, 1) - 127 + 7, 127);
    // output slots 4 lane .. 4 lane + 3 of the group, in MMA order
    uint32_t out[2] = {0, 0};
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        const int o = 4 * lane + j;
        int src, p;
        if (grid == kInt3) {
            const int ob = o & 31, r = ob >> 2, sl = ob & 3;
            const int f = kMmaFieldInt3[r][sl >> 1];
            src = (o & ~31) + 2 * f + (sl & 1);
            p = kPosInt3[f];
        } else {
            src = o;
            p = pos_int2((o & 15) >> 1);
        }
        const int sh = 133 - S - p;  // 1 .. 252: applied as two exact power-of-two factors
        const int s1 = sh >> 1, s2 = sh - s1;
        const float v = bf16_bits_to_float(xg[src]) * __int_as_float((s1 + 127) << 23) *
                        __int_as_float((s2 + 127) << 23);
        const uint32_t b = __bfloat16_as_ushort(__float2bfloat16_rn(v));  // exact: 8 significant bits
        out[j >> 1] |= b << (16 * (j & 1));
    }
    const float off = grid == kInt3 ? 4.f : 2.f;
    if (I.rec) {  // batch-1 record (M == 1)
        uint8_t* rec = I.rec + grp * kRecBytes;
        *reinterpret_cast<uint2*>(rec + 8 * lane + (lane >= 16 ? 16 : 0)) = make_uint2(out[0], out[1]);
        if (lane == 0)
            *reinterpret_cast<float4*>(rec + 128) = make_float4(off * sum, __int_as_float((S + 127) << 23), 0.f, 0.f);
        return;
    }
    *reinterpret_cast<uint2*>(I.xs + (int64_t)m * K + grp * kGroup + 4 * lane) = make_uint2(out[0], out[1]);
    if (lane == 0) I.cf[grp * M + m] = make_float2(off * sum, __int_as_float((S + 127) << 23));
}

// ---------------------------------------------------------------------------
// Main kernel.
//
// A warp owns a 32-row tile (two 16-row MMA tiles sharing every activation
// fragment) and a contiguous range of 128-groups of K; the item's ksplit (S)
// warps of a tile cover K and reduce in shared memory.  Shared memory per
// CTA: a ring of kStages group stages per warp (32 rows x one group of
// packed codes: 1 KB for 2 bits, 1.5 KB for 3), the warp's scales for its
// whole group range, and the cross-warp reduction buffer.
constexpr int kStages = 4;
constexpr int kStageBytes = 1536;
constexpr int kRingBytes = kWarps * kStages * kStageBytes;
constexpr int kRows = 32;  // rows per warp tile

template <int NT>
struct Cols {
    const uint16_t* xs[NT];   // prepared activations of column 8 nt + g, at 32 t of group gb
    const float2* cf[NT][2];  // (offset * sum, 2^S) of columns 8 nt + 2t, + 1, at group gb
};

template <int NT>
__device__ __forceinline__ void mma_tiles(float (&d)[2][NT][4], const uint32_t (&a)[2][4], const uint4 (&xv)[NT],
                                          bool hi) {
#pragma unroll
    for (int rt = 0; rt < 2; ++rt)
#pragma unroll
        for (int nt = 0; nt < NT; ++nt)
            mma16816(d[rt][nt], a[rt][0], a[rt][1], a[rt][2], a[rt][3], hi ? xv[nt].z : xv[nt].x,
                     hi ? xv[nt].w : xv[nt].y);
}

// One 128-group: decode the lane's codes of rows g, g+8 (MMA tile 0) and
// g+16, g+24 (MMA tile 1) from the stage, run the MMAs, scale, accumulate.
template <int KIND, int NT, bool M1>
__device__ __forceinline__ void group_step(const uint8_t* stage, int g, int t, const uint16_t* const (&xs)[NT],
                                           const float2* const (&cf)[NT][2], const float (&sc)[4],
                                           float (&acc)[2][NT][4]) {
    float d[2][NT][4];
#pragma unroll
    for (int rt = 0; rt < 2; ++rt)
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) d[rt][nt][0] = d[rt][nt][1] = d[rt][nt][2] = d[rt][nt][3] = 0.f;
    if (KIND == 0) {
        uint2 wv[4];
#pragma unroll
        for (int q = 0; q < 4; ++q) wv[q] = *reinterpret_cast<const uint2*>(stage + (g + 8 * q) * 32 + 8 * t);
#pragma unroll
        for (int w = 0; w < 2; ++w) {
            uint4 xv[2][NT];
#pragma unroll
            for (int nt = 0; nt < NT; ++nt) {
                xv[0][nt] = ld_act_u4(xs[nt] + 16 * w);
                xv[1][nt] = ld_act_u4(xs[nt] + 16 * w + 8);
            }
            uint32_t W[4], H[4];
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                W[q] = w ? wv[q].y : wv[q].x;
                H[q] = shr_fma(W[q], 8);
            }
#pragma unroll
            for (int r = 0; r < 4; ++r) {
                // fields 2r, 2r+1: r < 2 in place, r >= 2 from the >> 8 copy
                const uint32_t m0 = 0x00030003u << (4 * (r & 1)), m1 = 0x000C000Cu << (4 * (r & 1));
                uint32_t a[2][4];
#pragma unroll
                for (int rt = 0; rt < 2; ++rt) {
                    const uint32_t A = r < 2 ? W[2 * rt] : H[2 * rt], B = r < 2 ? W[2 * rt + 1] : H[2 * rt + 1];
                    a[rt][0] = A & m0;
                    a[rt][1] = B & m0;
                    a[rt][2] = A & m1;
                    a[rt][3] = B & m1;
                }
                mma_tiles<NT>(d, a, xv[r >> 1], r & 1);
            }
        }
    } else {
        uint32_t P[4][3];
#pragma unroll
        for (int q = 0; q < 4; ++q)
#pragma unroll
            for (int p = 0; p < 3; ++p)
                P[q][p] = *reinterpret_cast<const uint32_t*>(stage + (g + 8 * q) * 48 + 12 * t + 4 * p);
        uint4 xv[4][NT];
#pragma unroll
        for (int nt = 0; nt < NT; ++nt)
#pragma unroll
            for (int q = 0; q < 4; ++q) xv[q][nt] = ld_act_u4(xs[nt] + 8 * q);
        // planes 1 and 2 shifted left by 1 and 2: field m's three bits at m, m+1, m+2
        uint32_t q1[4], q2[4];
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            q1[q] = P[q][1] << 1;
            q2[q] = P[q][2] << 2;
        }
        uint32_t zA[4], zB[4];
#pragma unroll
        for (int q = 0; q < 4; ++q) {  // sets A (fields 0,3,6,9,12) and B (1,4,7,10,13)
            zA[q] = bit_mux(bit_mux(P[q][0], q1[q], bits_at(0, 5, 1)), q2[q], bits_at(0, 5, 2));
            zB[q] = bit_mux(bit_mux(P[q][0], q1[q], bits_at(1, 5, 1)), q2[q], bits_at(1, 5, 2));
        }
        auto emit = [&](int r, const uint32_t (&fa)[4], uint32_t ma, const uint32_t (&fb)[4], uint32_t mb) {
            uint32_t a[2][4];
#pragma unroll
            for (int rt = 0; rt < 2; ++rt) {
                a[rt][0] = fa[2 * rt] & ma;
                a[rt][1] = fa[2 * rt + 1] & ma;
                a[rt][2] = fb[2 * rt] & mb;
                a[rt][3] = fb[2 * rt + 1] & mb;
            }
            mma_tiles<NT>(d, a, xv[r >> 1], r & 1);
        };
        emit(0, zA, 0x00070007u, zB, 0x000E000Eu);
        emit(1, zA, 0x00380038u, zB, 0x00700070u);
        uint32_t s6A[4], s6B[4];
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            s6A[q] = shr_fma(zA[q], 6);
            s6B[q] = shr_fma(zB[q], 6);
        }
        emit(2, s6A, 0x00070007u, s6B, 0x000E000Eu);
        emit(3, s6A, 0x00380038u, s6B, 0x00700070u);
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            s6A[q] = shr_fma(zA[q], 12);
            s6B[q] = shr_fma(zB[q], 12);
        }
        emit(4, s6A, 0x00070007u, s6B, 0x000E000Eu);
        uint32_t zC[4], zC6[4];
#pragma unroll
        for (int q = 0; q < 4; ++q) {  // set C (fields 2,5,8,11)
            zC[q] = bit_mux(bit_mux(P[q][0], q1[q], bits_at(2, 4, 1)), q2[q], bits_at(2, 4, 2));
            zC6[q] = shr_fma(zC[q], 6);
        }
        emit(5, zC, 0x001C001Cu, zC, 0x00E000E0u);
        emit(6, zC6, 0x001C001Cu, zC6, 0x00E000E0u);
        // fields 14, 15 use plane bits 14/15 and 30/31, which the left shifts push out of the word:
        // realign the raw planes to the right instead, plane p by 14 - p, so plane p of field 14
        // lands at bit p (and 16 + p), of field 15 at bit p + 1 (and 17 + p)
        uint32_t z14[4], z15[4];
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            const uint32_t r0 = shr_fma(P[q][0], 14), r1 = shr_fma(P[q][1], 13), r2 = shr_fma(P[q][2], 12);
            z14[q] = bit_mux(bit_mux(r0, r1, 0x00020002u), r2, 0x00040004u);
            z15[q] = bit_mux(bit_mux(r0, r1, 0x00040004u), r2, 0x00080008u);
        }
        emit(7, z14, 0x00070007u, z15, 0x000E000Eu);
    }
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
        const float2 c0 = ld_act_f2(cf[nt][0]);
        const float2 c1 = M1 ? c0 : ld_act_f2(cf[nt][1]);
#pragma unroll
        for (int rt = 0; rt < 2; ++rt) {
            acc[rt][nt][0] = fmaf(sc[2 * rt], fmaf(c0.y, d[rt][nt][0], -c0.x), acc[rt][nt][0]);
            acc[rt][nt][2] = fmaf(sc[2 * rt + 1], fmaf(c0.y, d[rt][nt][2], -c0.x), acc[rt][nt][2]);
            if (!M1) {
                acc[rt][nt][1] = fmaf(sc[2 * rt], fmaf(c1.y, d[rt][nt][1], -c1.x), acc[rt][nt][1]);
                acc[rt][nt][3] = fmaf(sc[2 * rt + 1], fmaf(c1.y, d[rt][nt][3], -c1.x), acc[rt][nt][3]);
            }
        }
    }
}

template <int KIND, int NT, bool M1>
__device__ __forceinline__ void run_tile(const Item& I, int64_t cta_local, int scl_stride, uint8_t* smem) {
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int g = lane >> 2, t = lane & 3;
    const int S = I.ksplit;
    const int tl = warp / S, ks = warp - tl * S;
    const int64_t N = I.N, K = I.K, G = K / kGroup;
    const int M = I.M;
    const int64_t row0 = (cta_local * (kWarps / S) + tl) * kRows;
    const bool active = row0 < N;
    constexpr int RB = KIND == 0 ? 32 : 48;  // bytes of one row in one group
    const int64_t rbytes = KIND == 0 ? K / 4 : 3 * K / 8;
    const int64_t gb = G * ks / S, ge = G * (ks + 1) / S;
    const int ng = active ? (int)(ge - gb) : 0;

    uint8_t* ring = smem + warp * (kStages * kStageBytes);
    uint16_t* scl = reinterpret_cast<uint16_t*>(smem + kRingBytes) + warp * kRows * scl_stride;
    float* red = reinterpret_cast<float*>(smem + kRingBytes + kWarps * kRows * scl_stride * 2);

    // --- copies: the stage is kRows rows x RB bytes = (2 or 3) 16-byte chunks per lane;
    //     chunk c = lane + 32 i goes to row c / (RB/16), part c % (RB/16)
    constexpr int NCH = KIND == 0 ? 2 : 3;
    const uint8_t* src[NCH];
    uint32_t dst[NCH];
#pragma unroll
    for (int i = 0; i < NCH; ++i) {
        const int c = lane + 32 * i, r = c / (RB / 16), part = c % (RB / 16);
        const int64_t row = min(row0 + r, N - 1);
        src[i] = I.packed + row * rbytes + gb * RB + 16 * part;
        dst[i] = r * RB + 16 * part;
    }
    const uint32_t ring_s = smem_u32(ring);
    int issued = 0;
    auto issue = [&]() {  // copies of the warp's next group into stage issued % kStages
        if (issued < ng) {
            const uint32_t st = ring_s + (issued & (kStages - 1)) * kStageBytes;
#pragma unroll
            for (int i = 0; i < NCH; ++i) cp_async16(st + dst[i], src[i] + (int64_t)issued * RB);
        }
        ++issued;
        cp_commit();
    };
#pragma unroll
    for (int j = 0; j < kStages - 1; ++j) issue();

    // --- this warp's scales, all groups of its range: lane r stages row r (row r, group j at
    //     scl[r * stride + j]; stride = 2 mod 4 keeps the 32 rows in distinct banks)
    {
        const uint16_t* sp = I.scales + min(row0 + lane, N - 1) * G + gb;
        for (int j = 0; j < ng; ++j) scl[lane * scl_stride + j] = ld_stream_u16(sp + j);
    }

    const uint16_t* xs[NT];
    const float2* cf[NT][2];
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
        const int colB = nt * 8 + g, c0 = nt * 8 + 2 * t;
        xs[nt] = I.xs + (int64_t)(colB < M ? colB : M - 1) * K + 32 * t + gb * kGroup;
        cf[nt][0] = I.cf + (c0 < M ? c0 : M - 1) + gb * M;
        cf[nt][1] = I.cf + (c0 + 1 < M ? c0 + 1 : M - 1) + gb * M;
    }
    float acc[2][NT][4];
#pragma unroll
    for (int rt = 0; rt < 2; ++rt)
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) acc[rt][nt][0] = acc[rt][nt][1] = acc[rt][nt][2] = acc[rt][nt][3] = 0.f;

    pdl_wait();  // prepared activations are ready past this point
#pragma unroll 1
    for (int j = 0; j < ng; ++j) {
        cp_wait<kStages - 2>();
        __syncwarp();  // every lane's copies of this stage (and the scales) are visible
        const uint8_t* stage = ring + (j & (kStages - 1)) * kStageBytes;
        float sc[4];
#pragma unroll
        for (int q = 0; q < 4; ++q) sc[q] = bf16_bits_to_float(scl[(g + 8 * q) * scl_stride + j]);
        issue();  // refills the stage read in step j - 1 (every lane is past it)
        group_step<KIND, NT, M1>(stage, g, t, xs, cf, sc, acc);
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
            xs[nt] += kGroup;
            cf[nt][0] += M;
            cf[nt][1] += M;
        }
    }
    cp_wait<0>();

    constexpr int NV = 2 * NT * 4;  // accumulators per lane
    if (S > 1) {
#pragma unroll
        for (int rt = 0; rt < 2; ++rt)
#pragma unroll
            for (int nt = 0; nt < NT; ++nt)
#pragma unroll
                for (int i = 0; i < 4; ++i) red[(warp * NV + (rt * NT + nt) * 4 + i) * 32 + lane] = acc[rt][nt][i];
        __syncthreads();
        if (ks != 0 || !active) return;
#pragma unroll
        for (int rt = 0; rt < 2; ++rt)
#pragma unroll
            for (int nt = 0; nt < NT; ++nt)
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    float v = acc[rt][nt][i];
                    for (int s2 = 1; s2 < S; ++s2) v += red[((warp + s2) * NV + (rt * NT + nt) * 4 + i) * 32 + lane];
                    acc[rt][nt][i] = v;
                }
    } else if (!active) {
        return;
    }
#pragma unroll
    for (int rt = 0; rt < 2; ++rt)
#pragma unroll
        for (int nt = 0; nt < NT; ++nt)
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const int64_t row = row0 + 16 * rt + g + ((i >> 1) ? 8 : 0);
                const int col = nt * 8 + 2 * t + (i & 1);
                if (row < N && col < M && (!M1 || col == 0)) {
                    const float v = acc[rt][nt][i];
                    if (I.ydt == kF32) static_cast<float*>(I.Y)[(int64_t)col * I.ldy + row] = v;
                    else static_cast<__nv_bfloat16*>(I.Y)[(int64_t)col * I.ldy + row] = __float2bfloat16_rn(v);
                }
            }
}

template <int NT, bool M1>
__global__ void __launch_bounds__(kThreads, NT == 1 ? 3 : 2) k_linear(const __grid_constant__ Launch L) {
    extern __shared__ __align__(16) uint8_t smem[];
    // Every CTA of this grid is resident once all have passed this point, so
    // a dependent launch (the next overlapped call) cannot starve it.
    pdl_trigger();
    const int u = blockIdx.x;
    int ii = 0;
    for (int i = 1; i < L.n_items; ++i)
        if (u >= L.it[i].cta_begin) ii = i;
    const Item& I = L.it[ii];
    if (I.grid == kInt3) run_tile<1, NT, M1>(I, u - I.cta_begin, L.scl_stride, smem);
    else run_tile<0, NT, M1>(I, u - I.cta_begin, L.scl_stride, smem);
}

// ---------------------------------------------------------------------------
// Batch-1 kernel (k_gemv_tma): stream-K over TMA-staged chunks.
//
// Persistent warps, one contiguous equal-cost range of chunks each
// (tb_partition.h), across tile and item boundaries, so the copy ring never
// drains at a tile boundary.  A tile whose K the warp covers entirely is
// written directly; a tile shared by several warps is combined by the last
// of them to finish (per-tile arrival counter), which adds the partial sums
// in warp order, so the result does not depend on timing.
//
// Reading 32 rows x 32 bytes per warp with per-lane 16-byte copies leaves
// each load instruction touching 32 cache lines for 16 to 32 bytes apiece:
// on B200 that access pattern tops out near 4.5 TB/s however it is issued
// from the SM.  Here lane 0 of each warp instead issues one 2-D tensor copy
// per chunk -- 32 rows x 128 bytes (four 2-bit groups, 128-byte swizzled) or
// 32 rows x 96 bytes (two 3-bit groups) -- plus one bulk copy of the chunk's
// prepared activation records, into a two-stage ring; both complete on the
// stage's mbarrier.  Per group, the warp decodes its two 16-row MMA tiles
// with LOP3 masks and runs sixteen mma.sync m16n8k16 (bf16, fp32 accumulate).
constexpr int kTMStageB = 6144;                // weights box (<= 4 KB) + records (<= 4 x 272 B)
constexpr int kTMRec = 4096;                   // offset of the records in a stage
constexpr int kTMWarpB = 2 * kTMStageB;        // two stages per warp
constexpr int kTMSmem = kWarps * kTMWarpB + 1024;  // + alignment slack (swizzled boxes need 1 KB alignment)
constexpr long long kTMWaitCycles = 4000000000LL;  // about 2 s

__device__ unsigned int g_tm_timeouts = 0;  // bounded waits of k_gemv_tma that gave up

__device__ __forceinline__ void tm_bar_init(uint32_t bar) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;" ::"r"(bar) : "memory");
}
__device__ __forceinline__ void tm_expect(uint32_t bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes) : "memory");
}
// all lanes wait; true when the phase completed, false (counted) after about kTMWaitCycles
__device__ __forceinline__ bool tm_wait(uint32_t bar, uint32_t parity) {
    const long long t0 = clock64();
    for (;;) {
        uint32_t done;
        asm volatile(
            "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n selp.u32 %0, 1, 0, p;\n}"
            : "=r"(done)
            : "r"(bar), "r"(parity)
            : "memory");
        if (done) return true;
        if (clock64() - t0 > kTMWaitCycles) {
            atomicAdd(&g_tm_timeouts, 1u);
            return false;
        }
    }
}
// 2-D tiled tensor copy (no multicast): box at (x bytes, y rows) of map -> dst
__device__ __forceinline__ void tm_load_box(uint32_t dst, const CUtensorMap* map, int x, int y, uint32_t bar) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];" ::"r"(
            dst),
        "l"(map), "r"(x), "r"(y), "r"(bar)
        : "memory");
}
// 1-D bulk copy (no multicast)
__device__ __forceinline__ void tm_load_bulk(uint32_t dst, const void* src, uint32_t bytes, uint32_t bar) {
    asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(dst),
                 "l"(src), "r"(bytes), "r"(bar)
                 : "memory");
}

// One group gi of a chunk held in stage: 32 rows x 128 codes, two 16-row MMA
// tiles.  Weights: 2-bit rows are 128 bytes, 128-byte swizzled
// (16-byte unit u of row r at unit u ^ (r & 7)); 3-bit rows are 96 bytes.
template <int KIND>
__device__ __forceinline__ void tm_step(const uint8_t* stage, int gi, uint32_t srow, int g, int t, float (&acc)[4]) {
    float d[2][4];
    bool first = true;  // the first MMA of each chain starts from zero
    auto mma = [&](int rt, uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3, uint32_t b0, uint32_t b1) {
        if (first) mma16816_z(d[rt], a0, a1, a2, a3, b0, b1);
        else mma16816(d[rt], a0, a1, a2, a3, b0, b1);
    };
    const uint8_t* rec = stage + kTMRec + gi * kRecBytes;
    auto xfrag = [&](int q) {  // B fragment: codes 32 t + 8 q .. + 7 of the group
        const int c = 4 * t + q;
        return *reinterpret_cast<const uint4*>(rec + 16 * c + (c >= 8 ? 16 : 0));
    };
    if (KIND == 0) {
        uint2 wv[4];
        // row g + 8 q, bytes 32 gi + 8 t .. + 7: 16-byte unit 2 gi + t / 2, swizzled by (g + 8 q) & 7 = g
        const int off = (((2 * gi + (t >> 1)) ^ g) << 4) + 8 * (t & 1);
#pragma unroll
        for (int q = 0; q < 4; ++q) wv[q] = *reinterpret_cast<const uint2*>(stage + (g + 8 * q) * 128 + off);
#pragma unroll
        for (int w = 0; w < 2; ++w) {
            const uint4 xv0 = xfrag(2 * w), xv1 = xfrag(2 * w + 1);
            uint32_t W[4], H[4];
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                W[q] = w ? wv[q].y : wv[q].x;
                H[q] = shr_fma(W[q], 8);
            }
#pragma unroll
            for (int r = 0; r < 4; ++r) {
                const uint32_t m0 = 0x00030003u << (4 * (r & 1)), m1 = 0x000C000Cu << (4 * (r & 1));
                const uint4 v = (r >> 1) ? xv1 : xv0;
#pragma unroll
                for (int rt = 0; rt < 2; ++rt) {
                    const uint32_t A = r < 2 ? W[2 * rt] : H[2 * rt], B = r < 2 ? W[2 * rt + 1] : H[2 * rt + 1];
                    mma(rt, A & m0, B & m0, A & m1, B & m1, (r & 1) ? v.z : v.x, (r & 1) ? v.w : v.y);
                }
                first = false;
            }
        }
    } else {
        uint4 xv[4];
#pragma unroll
        for (int q = 0; q < 4; ++q) xv[q] = xfrag(q);
#pragma unroll
        for (int rt = 0; rt < 2; ++rt) {
            uint32_t P[2][3];
#pragma unroll
            for (int h = 0; h < 2; ++h)
#pragma unroll
                for (int p = 0; p < 3; ++p)
                    P[h][p] = *reinterpret_cast<const uint32_t*>(stage + (g + 8 * (2 * rt + h)) * 96 + 48 * gi + 12 * t +
                                                                 4 * p);
            uint32_t q1[2], q2[2], zA[2], zB[2];
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                q1[h] = P[h][1] << 1;
                q2[h] = P[h][2] << 2;
                zA[h] = bit_mux(bit_mux(P[h][0], q1[h], bits_at(0, 5, 1)), q2[h], bits_at(0, 5, 2));
                zB[h] = bit_mux(bit_mux(P[h][0], q1[h], bits_at(1, 5, 1)), q2[h], bits_at(1, 5, 2));
            }
            bool first3 = true;
            auto emit = [&](int r, const uint32_t (&fa)[2], uint32_t ma, const uint32_t (&fb)[2], uint32_t mb) {
                const uint4 v = xv[r >> 1];
                if (first3) mma16816_z(d[rt], fa[0] & ma, fa[1] & ma, fb[0] & mb, fb[1] & mb, (r & 1) ? v.z : v.x,
                                       (r & 1) ? v.w : v.y);
                else mma16816(d[rt], fa[0] & ma, fa[1] & ma, fb[0] & mb, fb[1] & mb, (r & 1) ? v.z : v.x,
                              (r & 1) ? v.w : v.y);
                first3 = false;
            };
            emit(0, zA, 0x00070007u, zB, 0x000E000Eu);
            emit(1, zA, 0x00380038u, zB, 0x00700070u);
            uint32_t sA[2], sB[2];
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                sA[h] = shr_fma(zA[h], 6);
                sB[h] = shr_fma(zB[h], 6);
            }
            emit(2, sA, 0x00070007u, sB, 0x000E000Eu);
            emit(3, sA, 0x00380038u, sB, 0x00700070u);
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                sA[h] = shr_fma(zA[h], 12);
                sB[h] = shr_fma(zB[h], 12);
            }
            emit(4, sA, 0x00070007u, sB, 0x000E000Eu);
            uint32_t zC[2], zC6[2];
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                zC[h] = bit_mux(bit_mux(P[h][0], q1[h], bits_at(2, 4, 1)), q2[h], bits_at(2, 4, 2));
                zC6[h] = shr_fma(zC[h], 6);
            }
            emit(5, zC, 0x001C001Cu, zC, 0x00E000E0u);
            emit(6, zC6, 0x001C001Cu, zC6, 0x00E000E0u);
            uint32_t z14[2], z15[2];
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                const uint32_t r0 = shr_fma(P[h][0], 14), r1 = shr_fma(P[h][1], 13), r2 = shr_fma(P[h][2], 12);
                z14[h] = bit_mux(bit_mux(r0, r1, 0x00020002u), r2, 0x00040004u);
                z15[h] = bit_mux(bit_mux(r0, r1, 0x00040004u), r2, 0x00080008u);
            }
            emit(7, z14, 0x00070007u, z15, 0x000E000Eu);
        }
    }
    const float2 c = *reinterpret_cast<const float2*>(rec + 128);
    float sc[4];
#pragma unroll
    for (int q = 0; q < 4; ++q) sc[q] = bf16_bits_to_float(__shfl_sync(0xffffffffu, srow, g + 8 * q));
#pragma unroll
    for (int rt = 0; rt < 2; ++rt) {
        acc[2 * rt] = fmaf(sc[2 * rt], fmaf(c.y, d[rt][0], -c.x), acc[2 * rt]);
        acc[2 * rt + 1] = fmaf(sc[2 * rt + 1], fmaf(c.y, d[rt][2], -c.x), acc[2 * rt + 1]);
    }
}

// End of a warp's segment of a tile: write y, or hand the partial sums over
// and combine them if this warp arrives last (the contributors
// are the owners of the tile's first and last chunk start -- every warp in
// between owns at least one chunk start because the launcher keeps the
// quota at least one chunk's cost).
__device__ __noinline__ void tm_flush(const TMLaunch& L, int part, int64_t wg, int item, uint32_t tile, bool whole,
                                      bool first_seg, float v0, float v1, float v2, float v3) {
    const TMItem& I = L.it[item];
    const SKPart& P = L.part[part];
    const int lane = threadIdx.x & 31, g = lane >> 2, t = lane & 3;
    const int64_t row0 = (int64_t)tile * kRows;
    const float v[4] = {v0, v1, v2, v3};
    if (whole) {
        if (t == 0) {
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                const int64_t row = row0 + g + 8 * q;
                if (row < I.N) {
                    if (I.ydt == kF32) static_cast<float*>(I.Y)[row] = v[q];
                    else static_cast<__nv_bfloat16*>(I.Y)[row] = __float2bfloat16_rn(v[q]);
                }
            }
        }
        return;
    }
    float* mine = L.partials + (wg * 2 + (first_seg ? 0 : 1)) * kRows;
    if (t == 0) {
#pragma unroll
        for (int q = 0; q < 4; ++q) __stcg(mine + g + 8 * q, v[q]);
    }
    __threadfence();
    __syncwarp();
    const uint32_t uc = (uint32_t)I.unit_cost;
    const uint32_t pA = (uint32_t)I.cost_base + tile * (uint32_t)I.G * uc;
    const uint32_t pZ = pA + (uint32_t)(I.cpt - 1) * (uint32_t)I.C * uc;
    const uint32_t w0 = part_owner(pA, P.Q), w1 = part_owner(pZ, P.Q);
    int last = 0;
    if (lane == 0) last = atomicAdd(L.counters + I.tile_base + tile, 1) == (int)(w1 - w0);
    last = __shfl_sync(0xffffffffu, last, 0);
    if (!last) return;
    __threadfence();
    const uint32_t cA = (uint32_t)I.chunk_base + tile * (uint32_t)I.cpt;
    float sum = 0.f;
    for (uint32_t w = w0; w <= w1; ++w) {
        // a warp that starts inside this tile has it as its first segment (slot 0), an earlier one
        // as its last (slot 1)
        const uint32_t wb = part_first_chunk(L.it + P.first, P.count, w * P.Q);
        sum += __ldcg(L.partials + ((int64_t)(P.W0 + w) * 2 + (wb >= cA ? 0 : 1)) * kRows + lane);
    }
    const int64_t row = row0 + lane;
    if (row < I.N) {
        if (I.ydt == kF32) static_cast<float*>(I.Y)[row] = sum;
        else static_cast<__nv_bfloat16*>(I.Y)[row] = __float2bfloat16_rn(sum);
    }
}

// One warp of k_gemv_tma for code width KIND (0: 2-bit container, 1: 3-bit).
template <int KIND>
__device__ __forceinline__ void tm_warp(const TMLaunch& L, int part, uint32_t w, int64_t wg, uint8_t* base,
                                        uint64_t* bars) {
    constexpr int C = KIND ? 2 : 4;         // groups per chunk
    constexpr int WB = C * (KIND ? 48 : 32);  // box width in bytes: 96 or 128
    const SKPart& P = L.part[part];
    const TMItem* items = L.it + P.first;
    const CUtensorMap* maps = L.maps + P.first;
    const int lane = threadIdx.x & 31, g = lane >> 2, t = lane & 3;
    uint32_t cb, ce;
    part_chunk_range(items, P.count, w, P.Q, P.C, &cb, &ce);
    if (cb >= ce) return;
    const int32_t n = (int32_t)(ce - cb);
    const uint32_t base_s = smem_u32(base);
    const uint32_t bar0 = smem_u32(bars), bar1 = bar0 + 8;

    // ---- locate the first chunk
    int c_item = 0;
    for (int i = 1; i < P.count; ++i)
        if (cb >= (uint32_t)items[i].chunk_base) c_item = i;
    uint32_t c_tile;
    int32_t c_j;
    {
        const uint32_t local = cb - (uint32_t)items[c_item].chunk_base, cpt = (uint32_t)items[c_item].cpt;
        c_tile = local / cpt;
        c_j = (int32_t)(local - c_tile * cpt);
    }

    // The fields of the item under each cursor live in registers and are
    // re-read (from the kernel parameters, through a dynamic index) only when
    // the cursor moves on to another item.
    struct Cur {
        const uint16_t* scales;
        const uint8_t* rec;
        int64_t N;
        int32_t G, cpt, T;
    };
    auto cur_of = [&](int i) {
        const TMItem& I = items[i];
        return Cur{I.scales, I.rec, I.N, I.G, I.cpt, I.T};
    };

    // ---- issue cursor: lane 0 copies, every lane loads its row's scales
    int i_item = c_item;
    uint32_t i_tile = c_tile;
    int32_t i_j = c_j;
    Cur ic = cur_of(i_item);
    auto issue = [&](uint32_t st, uint32_t bar, bool box, bool recs, uint32_t (&sc)[C]) {
        const int geff = min(C, ic.G - i_j * C);
        if (lane == 0) {
            if (box) {
                asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
                tm_expect(bar, (uint32_t)(32 * WB + geff * kRecBytes));
                tm_load_box(st, &maps[i_item], i_j * WB, (int)(i_tile * kRows), bar);
            }
            if (recs) tm_load_bulk(st + kTMRec, ic.rec + (int64_t)i_j * C * kRecBytes, (uint32_t)(geff * kRecBytes), bar);
        }
        if (box) {
            const int64_t row = min((int64_t)i_tile * kRows + lane, ic.N - 1);
            const uint16_t* sp = ic.scales + row * ic.G + i_j * C;
#pragma unroll
            for (int k = 0; k < C; ++k) sc[k] = k < geff ? (uint32_t)__ldg(sp + k) : 0u;
        }
    };
    auto advance = [&]() {
        if (++i_j == ic.cpt) {
            i_j = 0;
            if (++i_tile == (uint32_t)ic.T) {
                i_tile = 0;
                if (++i_item < P.count) ic = cur_of(i_item);
            }
        }
    };

    uint32_t sc[2][C];
    // first chunk: weights and scales before the preparation kernel is waited for, records after
    issue(base_s, bar0, true, false, sc[0]);
    pdl_wait();  // prepared records and zeroed tile counters are ready past this point
    issue(base_s, bar0, false, true, sc[0]);
    advance();

    int32_t seg_j = c_j;
    bool first_seg = true;
    Cur cc = cur_of(c_item);
    float acc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll 1
    for (int32_t k0 = 0; k0 < n; k0 += 2) {
#pragma unroll
        for (int u = 0; u < 2; ++u) {
            const int32_t k = k0 + u;
            if (k < n) {
                // stage 1 - u held chunk k - 1, which every lane finished (syncwarp below)
                if (k + 1 < n) {
                    issue(base_s + (1 - u) * kTMStageB, u ? bar0 : bar1, true, true, sc[1 - u]);
                    advance();
                }
                if (!__all_sync(0xffffffffu, tm_wait(u ? bar1 : bar0, (uint32_t)(k >> 1) & 1u))) {
                    // give up: let the other stage's copy land (bounded) before leaving
                    if (k + 1 < n) tm_wait(u ? bar0 : bar1, (uint32_t)((k + 1) >> 1) & 1u);
                    return;
                }
                const uint8_t* stage = base + u * kTMStageB;
                const int geff = min(C, cc.G - c_j * C);
#pragma unroll
                for (int gi = 0; gi < C; ++gi)
                    if (gi < geff) tm_step<KIND>(stage, gi, sc[u][gi], g, t, acc);
                ++c_j;
                const bool more = k + 1 < n;
                if (c_j == cc.cpt || !more) {
                    tm_flush(L, part, wg, P.first + c_item, c_tile, seg_j == 0 && c_j == cc.cpt, first_seg, acc[0],
                             acc[1], acc[2], acc[3]);
                    acc[0] = acc[1] = acc[2] = acc[3] = 0.f;
                    first_seg = false;
                    seg_j = c_j = 0;
                    if (more && ++c_tile == (uint32_t)cc.T) {
                        c_tile = 0;
                        cc = cur_of(++c_item);  // more chunks follow, so the next item exists
                    }
                }
                __syncwarp();
            }
        }
    }
}

__global__ void __launch_bounds__(kThreads, 2) k_gemv_tma(const __grid_constant__ TMLaunch L) {
    extern __shared__ uint8_t smem_raw[];
    __shared__ __align__(8) uint64_t bars[kWarps][2];
    pdl_trigger();
    const int warp = threadIdx.x >> 5;
    const int64_t wg = (int64_t)blockIdx.x * kWarps + warp;
    if (wg >= L.W) return;  // whole warps; the kernel has no CTA-wide barrier
    // stages start on 1 KB boundaries (the 128-byte swizzle pattern repeats every 1 KB)
    const uint32_t raw = smem_u32(smem_raw);
    uint8_t* base = smem_raw + (((raw + 1023u) & ~1023u) - raw) + warp * kTMWarpB;
    if ((threadIdx.x & 31) == 0) {
        tm_bar_init(smem_u32(&bars[warp][0]));
        tm_bar_init(smem_u32(&bars[warp][1]));
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    __syncwarp();
    if (wg < L.part[0].W0 + L.part[0].W) tm_warp<1>(L, 0, (uint32_t)(wg - L.part[0].W0), wg, base, bars[warp]);
    else tm_warp<0>(L, 1, (uint32_t)(wg - L.part[1].W0), wg, base, bars[warp]);
}

cudaError_t launch_pdl(const void* fn, void** args, unsigned grid, size_t smem, cudaStream_t st, bool pdl) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(grid);
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = pdl ? 1 : 0;
    return cudaLaunchKernelExC(&cfg, fn, args);
}

// The dynamic shared memory limit is raised once per device and kernel (to
// the largest size any launch may ask for), so that later launches, including
// ones recorded into a CUDA graph, make no attribute calls.
template <int NT, bool M1>
cudaError_t launch_main(const Launch& L, int ctas, size_t smem, cudaStream_t st) {
    const void* fn = (const void*)k_linear<NT, M1>;
    static bool ready[64] = {false};
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= 64 || !ready[dev]) {
        e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, 227 * 1024);
        if (e != cudaSuccess) return e;
        if (dev >= 0 && dev < 64) ready[dev] = true;
    }
    void* args[] = {const_cast<Launch*>(&L)};
    return launch_pdl(fn, args, (unsigned)ctas, smem, st, true);
}


// ---- batch-1 TMA kernel: host side -------------------------------------------

typedef CUresult (*TMEncodeFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                               const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                               CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

// the driver's tensor-map encoder, looked up once through the runtime
TMEncodeFn tm_encoder() {
    static TMEncodeFn fn = []() -> TMEncodeFn {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) != cudaSuccess ||
            q != cudaDriverEntryPointSuccess)
            return nullptr;
        return reinterpret_cast<TMEncodeFn>(p);
    }();
    return fn;
}

bool tm_prepare_device(int dev) {
    static bool ready[64] = {false};
    if (dev < 0 || dev >= 64) return false;
    if (!ready[dev]) {
        if (cudaFuncSetAttribute((const void*)k_gemv_tma, cudaFuncAttributeMaxDynamicSharedMemorySize, kTMSmem) !=
            cudaSuccess)
            return false;
        ready[dev] = true;
    }
    return true;
}

}  // namespace

// Tensor map of one packed matrix for k_gemv_tma: bytes x rows, box of one
// chunk (128 bytes = four 2-bit groups, 128-byte swizzled; 96 bytes = two
// 3-bit groups) x 32 rows; rows and bytes past the end read as zero.
bool encode_gemv_tma_map(CUtensorMap* map, const void* packed, int grid, int64_t N, int64_t K) {
    TMEncodeFn enc = tm_encoder();
    if (!enc) return false;
    const bool three = grid == kInt3;
    const cuuint64_t dims[2] = {(cuuint64_t)row_bytes(grid, K), (cuuint64_t)N};
    const cuuint64_t strides[1] = {(cuuint64_t)row_bytes(grid, K)};
    const cuuint32_t box[2] = {three ? 96u : 128u, (cuuint32_t)kRows};
    const cuuint32_t es[2] = {1, 1};
    return enc(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(packed), dims, strides, box, es,
               CU_TENSOR_MAP_INTERLEAVE_NONE, three ? CU_TENSOR_MAP_SWIZZLE_NONE : CU_TENSOR_MAP_SWIZZLE_128B,
               CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

cudaError_t launch_gemv_tma(const Launch& P, int prep_warps, const TMLaunch& L, int ctas, bool overlap,
                            cudaStream_t st) {
    {
        void* args[] = {const_cast<Launch*>(&P), &prep_warps};
        cudaError_t e = launch_pdl((const void*)k_prep, args,
                                   (unsigned)std::max((prep_warps + kWarps - 1) / kWarps, 1), 0, st, overlap);
        if (e != cudaSuccess) return e;
    }
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (!tm_prepare_device(dev)) return cudaErrorInvalidDevice;
    void* args[] = {const_cast<TMLaunch*>(&L)};
    return launch_pdl((const void*)k_gemv_tma, args, (unsigned)ctas, kTMSmem, st, true);
}

// Warps of k_gemv_tma resident at once on the current device.
int gemv_tma_resident_warps() {
    static int warps[64] = {0};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 0;
    if (warps[dev] == 0) {
        int sms = 0, per_sm = 0;
        if (!tm_prepare_device(dev)) return 0;
        if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return 0;
        if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, k_gemv_tma, kThreads, kTMSmem) != cudaSuccess ||
            per_sm < 1)
            return 0;
        warps[dev] = sms * per_sm * kWarps;
    }
    return warps[dev];
}

unsigned int take_gemv_timeouts() {
    unsigned int v = 0, z = 0;
    if (cudaMemcpyFromSymbol(&v, g_tm_timeouts, sizeof(v)) != cudaSuccess) return 0xFFFFFFFFu;
    if (cudaMemcpyToSymbol(g_tm_timeouts, &z, sizeof(z)) != cudaSuccess) return 0xFFFFFFFFu;
    return v;
}

size_t linear_smem_bytes(int nt, int scl_stride) {
    return (size_t)kRingBytes + (size_t)kWarps * kRows * scl_stride * 2 + (size_t)kWarps * 2 * nt * 4 * 32 * 4;
}

cudaError_t launch_linear(const Launch& L, int nt, int ctas, int prep_warps, bool overlap, cudaStream_t st) {
    {
        void* args[] = {const_cast<Launch*>(&L), &prep_warps};
        cudaError_t e = launch_pdl((const void*)k_prep, args, (unsigned)((prep_warps + kWarps - 1) / kWarps), 0,
                                   st, overlap);
        if (e != cudaSuccess) return e;
    }
    bool m1 = true;
    for (int i = 0; i < L.n_items; ++i) m1 = m1 && L.it[i].M == 1;
    const size_t smem = linear_smem_bytes(nt, L.scl_stride);
    if (nt == 1) return m1 ? launch_main<1, true>(L, ctas, smem, st) : launch_main<1, false>(L, ctas, smem, st);
    return launch_main<2, false>(L, ctas, smem, st);
}

}  // namespace tb
