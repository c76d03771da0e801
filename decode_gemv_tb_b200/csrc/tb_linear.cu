// tb_linear.cu -- Y = X W^T for small batches (2 <= M <= 16 rows per
// launch) straight from the packed 2- and 3-bit codewords.
//
// ThinkBit page "ThinkBit은 2비트 양자화에서 추론 능력 보존을 추론 평가로
// 검증한다" (onedev.kr/papers/1416): section 어떻게 동작하나 -- w = c * s, one
// bf16 scale per 128 weights, dequantization is one multiply; section
// 무엇인가 -- decode reads every weight, so at small batch the product is
// bound by memory bandwidth.
//
// The arithmetic per output row n, batch row m and 128-group g is
//     Y[m][n] += s[n][g] * sum_k c[n][k] X[m][k]
// with the codeword c decoded exactly to bf16 (tb_device.cuh: the stored
// field OR'ed into the mantissa of 2^(7-p), minus 2^(7-p) + offset, two
// codes per LOP3 and one bf16x2 subtraction), so the tensor cores (mma.sync
// m16n8k16, bf16 in, fp32 accumulate) form every product c * x exactly and a
// zero codeword contributes nothing.  The decode keeps the codes in their
// natural order, so the B fragments are the activations themselves, read
// from X as they are (no preparation kernel, no workspace).
//
// Work split: a CTA of 8 warps owns 8/S tiles of 32 rows; the S warps of a
// tile split K by contiguous 128-groups and reduce through shared memory in
// a fixed order (deterministic, no atomics).  Each warp streams its rows'
// packed codes into a private shared-memory ring with L1-bypassing cp.async
// copies, kStages - 1 groups ahead.
#include "tb_device.cuh"
#include "tb_internal.h"

#include <algorithm>

namespace tb {
namespace {

constexpr int kWarps = 8;
constexpr int kThreads = kWarps * 32;

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
// A warp owns a 32-row tile (two 16-row MMA tiles sharing every activation
// fragment) and a contiguous range of 128-groups of K; the item's ksplit (S)
// warps of a tile cover K and reduce in shared memory.  Shared memory per
// CTA: a ring of kStages group stages per warp (32 rows x one group of
// packed codes: 1 KB for 2 bits, 1.5 KB for 3), the warp's scales for its
// whole group range, and the cross-warp reduction buffer.
//
// Lane (g, t) decodes codes 32t .. 32t+31 of each group of rows g, g+8
// (MMA tile 0) and g+16, g+24 (tile 1): two 2-bit words or one 3-bit plane
// triple per row, as sixteen bf16 pairs in natural order.  MMA i (0..7)
// takes pair 2i (codes 32t+4i, +1) in k slots 2t, 2t+1 and pair 2i+1
// (codes 32t+4i+2, +3) in slots 2t+8, 2t+9, so its B fragment is
// X[m][32t+4i .. 32t+4i+3]: the lane reads X[m][32t .. 32t+31] of the group,
// 64 contiguous bytes.
constexpr int kStages = 4;
constexpr int kStageBytes = 1536;
constexpr int kRingBytes = kWarps * kStages * kStageBytes;
constexpr int kRows = 32;  // rows per warp tile

template <int NT>
__device__ __forceinline__ void mma_pairs(float (&d)[2][NT][4], const uint32_t (&a)[2][4], const uint4 (&xv)[NT],
                                          bool hi) {
#pragma unroll
    for (int rt = 0; rt < 2; ++rt)
#pragma unroll
        for (int nt = 0; nt < NT; ++nt)
            mma16816(d[rt][nt], a[rt][0], a[rt][1], a[rt][2], a[rt][3], hi ? xv[nt].z : xv[nt].x,
                     hi ? xv[nt].w : xv[nt].y);
}

// One 128-group: decode the lane's codes of its four rows from the stage,
// run the MMAs, scale, accumulate.
template <int KIND, int NT>
__device__ __forceinline__ void group_step(const uint8_t* stage, int g, int t, const uint16_t* const (&xg)[NT],
                                           const float (&sc)[4], float (&acc)[2][NT][4]) {
    float d[2][NT][4];
#pragma unroll
    for (int rt = 0; rt < 2; ++rt)
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) d[rt][nt][0] = d[rt][nt][1] = d[rt][nt][2] = d[rt][nt][3] = 0.f;
    if (KIND == 0) {
        uint2 wv[4];  // row g + 8 q: words 2t, 2t+1 of the group
#pragma unroll
        for (int q = 0; q < 4; ++q) wv[q] = *reinterpret_cast<const uint2*>(stage + (g + 8 * q) * 32 + 8 * t);
#pragma unroll
        for (int w = 0; w < 2; ++w) {  // word w: codes 32t + 16w .. + 15, MMAs 4w .. 4w+3
            uint32_t r[4][8];
#pragma unroll
            for (int q = 0; q < 4; ++q) decode2_signed<2>(w ? wv[q].y : wv[q].x, r[q]);
#pragma unroll
            for (int h = 0; h < 2; ++h) {  // x[32t + 16w + 8h .. + 7]: MMAs 4w + 2h, 4w + 2h + 1
                uint4 xv[NT];
#pragma unroll
                for (int nt = 0; nt < NT; ++nt) xv[nt] = ld_act_u4(xg[nt] + 16 * w + 8 * h);
#pragma unroll
                for (int e = 0; e < 2; ++e) {
                    const int f = 4 * h + 2 * e;  // pairs f, f+1 of the word
                    const uint32_t a[2][4] = {{r[0][f], r[1][f], r[0][f + 1], r[1][f + 1]},
                                              {r[2][f], r[3][f], r[2][f + 1], r[3][f + 1]}};
                    mma_pairs<NT>(d, a, xv, e != 0);
                }
            }
        }
    } else {
        uint32_t r[4][16];  // row g + 8 q: the plane triple at bytes 12t of the group
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            const uint32_t* p = reinterpret_cast<const uint32_t*>(stage + (g + 8 * q) * 48 + 12 * t);
            decode3_signed(p[0], p[1], p[2], r[q]);
        }
#pragma unroll
        for (int h = 0; h < 4; ++h) {  // x[32t + 8h .. + 7]: MMAs 2h, 2h + 1
            uint4 xv[NT];
#pragma unroll
            for (int nt = 0; nt < NT; ++nt) xv[nt] = ld_act_u4(xg[nt] + 8 * h);
#pragma unroll
            for (int e = 0; e < 2; ++e) {
                const int f = 4 * h + 2 * e;
                const uint32_t a[2][4] = {{r[0][f], r[1][f], r[0][f + 1], r[1][f + 1]},
                                          {r[2][f], r[3][f], r[2][f + 1], r[3][f + 1]}};
                mma_pairs<NT>(d, a, xv, e != 0);
            }
        }
    }
#pragma unroll
    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
        for (int rt = 0; rt < 2; ++rt) {
            acc[rt][nt][0] = fmaf(sc[2 * rt], d[rt][nt][0], acc[rt][nt][0]);
            acc[rt][nt][1] = fmaf(sc[2 * rt], d[rt][nt][1], acc[rt][nt][1]);
            acc[rt][nt][2] = fmaf(sc[2 * rt + 1], d[rt][nt][2], acc[rt][nt][2]);
            acc[rt][nt][3] = fmaf(sc[2 * rt + 1], d[rt][nt][3], acc[rt][nt][3]);
        }
}

template <int KIND, int NT>
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

    // activations of batch row 8 nt + g (clamped: rows past M are computed and dropped)
    const uint16_t* xg[NT];
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
        const int m = nt * 8 + g;
        xg[nt] = I.X + (int64_t)(m < M ? m : M - 1) * I.ldx + gb * kGroup + 32 * t;
    }
    float acc[2][NT][4];
#pragma unroll
    for (int rt = 0; rt < 2; ++rt)
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) acc[rt][nt][0] = acc[rt][nt][1] = acc[rt][nt][2] = acc[rt][nt][3] = 0.f;

#pragma unroll 1
    for (int j = 0; j < ng; ++j) {
        cp_wait<kStages - 2>();
        __syncwarp();  // every lane's copies of this stage (and the scales) are visible
        const uint8_t* stage = ring + (j & (kStages - 1)) * kStageBytes;
        float sc[4];
#pragma unroll
        for (int q = 0; q < 4; ++q) sc[q] = bf16_bits_to_float(scl[(g + 8 * q) * scl_stride + j]);
        issue();  // refills the stage read in step j - 1 (every lane is past it)
        group_step<KIND, NT>(stage, g, t, xg, sc, acc);
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) xg[nt] += kGroup;
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
                if (row < N && col < M) {
                    const float v = acc[rt][nt][i];
                    if (I.ydt == kF32) static_cast<float*>(I.Y)[(int64_t)col * I.ldy + row] = v;
                    else static_cast<__nv_bfloat16*>(I.Y)[(int64_t)col * I.ldy + row] = __float2bfloat16_rn(v);
                }
            }
}

template <int NT>
__global__ void __launch_bounds__(kThreads, 2) k_linear(const __grid_constant__ Launch L) {
    extern __shared__ __align__(16) uint8_t smem[];
    const int u = blockIdx.x;
    int ii = 0;
    for (int i = 1; i < L.n_items; ++i)
        if (u >= L.it[i].cta_begin) ii = i;
    const Item& I = L.it[ii];
    if (I.grid == kInt3) run_tile<1, NT>(I, u - I.cta_begin, L.scl_stride, smem);
    else run_tile<0, NT>(I, u - I.cta_begin, L.scl_stride, smem);
}

// The dynamic shared memory limit is raised once per device and kernel (to
// the largest size any launch may ask for), so that later launches, including
// ones recorded into a CUDA graph, make no attribute calls.
template <int NT>
cudaError_t launch_main(const Launch& L, int ctas, size_t smem, cudaStream_t st) {
    const void* fn = (const void*)k_linear<NT>;
    static bool ready[64] = {false};
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= 64 || !ready[dev]) {
        e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, 227 * 1024);
        if (e != cudaSuccess) return e;
        if (dev >= 0 && dev < 64) ready[dev] = true;
    }
    k_linear<NT><<<(unsigned)ctas, kThreads, smem, st>>>(L);
    return cudaGetLastError();
}

}  // namespace

size_t linear_smem_bytes(int nt, int scl_stride) {
    return (size_t)kRingBytes + (size_t)kWarps * kRows * scl_stride * 2 + (size_t)kWarps * 2 * nt * 4 * 32 * 4;
}

cudaError_t launch_linear(const Launch& L, int nt, int ctas, cudaStream_t st) {
    const size_t smem = linear_smem_bytes(nt, L.scl_stride);
    return nt == 1 ? launch_main<1>(L, ctas, smem, st) : launch_main<2>(L, ctas, smem, st);
}

}  // namespace tb
