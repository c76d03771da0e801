// tb_pack.cu -- group scales, round-to-nearest quantize + bit-pack, unpack.
//
// ThinkBit page "ThinkBit은 2비트 양자화에서 추론 능력 보존을 추론 평가로
// 검증한다" (onedev.kr/papers/1416), section 어떻게 동작하나: w = c * s with
// one bf16 scale per 128 weights and a per-layer grid; section 무엇과
// 다른가: codewords are produced by rounding.  Tie rule, scale rule and the
// bit layout are the library's (include/tb.h).
//
// The 5-trits-per-byte ternary layout has its own pack and unpack kernels.
// All of them are HBM-bound streams: scales read the weights once,
// pack reads weights + scales and writes the packed codes, unpack reads
// the codes and writes one int8 per weight.
#include "tb_device.cuh"
#include "tb_internal.h"

namespace tb {
namespace {

// ---- weight loads -----------------------------------------------------------
template <int WT>
struct WLoad;
template <>
struct WLoad<kF32> {
    // 4 consecutive fp32
    static __device__ __forceinline__ void four(const void* base, int64_t idx, float (&v)[4]) {
        float4 f = __ldg(reinterpret_cast<const float4*>(static_cast<const float*>(base) + idx));
        v[0] = f.x; v[1] = f.y; v[2] = f.z; v[3] = f.w;
    }
    static __device__ __forceinline__ float one(const void* base, int64_t idx) {
        return __ldg(static_cast<const float*>(base) + idx);
    }
};
template <>
struct WLoad<kBF16> {
    static __device__ __forceinline__ void four(const void* base, int64_t idx, float (&v)[4]) {
        uint2 h = __ldg(reinterpret_cast<const uint2*>(static_cast<const uint16_t*>(base) + idx));
        v[0] = __uint_as_float(h.x << 16);
        v[1] = __uint_as_float(h.x & 0xFFFF0000u);
        v[2] = __uint_as_float(h.y << 16);
        v[3] = __uint_as_float(h.y & 0xFFFF0000u);
    }
    static __device__ __forceinline__ float one(const void* base, int64_t idx) {
        return __uint_as_float((uint32_t)__ldg(static_cast<const uint16_t*>(base) + idx) << 16);
    }
};

// ---- scales: one warp per (row, group) ---------------------------------------
template <int WT>
__global__ void __launch_bounds__(256) k_scales(const void* __restrict__ W, int64_t N, int64_t K, int grid,
                                                uint16_t* __restrict__ S) {
    const int64_t G = K / kGroup;
    const int64_t gw = (int64_t)blockIdx.x * 8 + (threadIdx.x >> 5);
    const int lane = threadIdx.x & 31;
    if (gw >= N * G) return;
    const int64_t n = gw / G, j = gw - n * G;
    float v[4];
    WLoad<WT>::four(W, n * K + j * kGroup + 4 * lane, v);
    float m = 0.f;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        float a = fabsf(v[i]);
        m = (a <= 3.402823466e38f) ? fmaxf(m, a) : m;  // finite entries only (NaN fails the compare)
    }
#pragma unroll
    for (int o = 16; o; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
    if (lane == 0) {
        // absmax / |qmin|, |qmin| a power of two: the product is the exact quotient, rounded once
        const float inv_d = grid == kTernary ? 1.f : (grid == kInt2 ? 0.5f : 0.25f);
        uint16_t s = __bfloat16_as_ushort(__float2bfloat16_rn(m * inv_d));
        if ((s & 0x7FFFu) == 0) s = 0x3F80;       // zero scale -> 1.0
        if ((s & 0x7FFFu) == 0x7F80u) s = 0x7F7F; // infinite scale -> largest finite bf16
        S[gw] = s;
    }
}

// ---- exact round-half-even quantization ------------------------------------------
// Per-group scale state.  mode 0: invalid scale (code 0, counted);
// mode 1: normal; mode 2: tiny scale, both operands pre-scaled by 2^64 so
// the residuals below never underflow.
struct QScale {
    float s, r;
    int mode;
};

__device__ __forceinline__ QScale make_qscale(uint16_t sbits) {
    QScale q;
    float s = bf16_bits_to_float(sbits);
    if (!(s > 0.f) || !(s <= 3.402823466e38f)) {
        q.mode = 0; q.s = 1.f; q.r = 1.f;
    } else if (s < 0x1p-60f) {
        q.mode = 2; q.s = s * 0x1p64f; q.r = 1.f / q.s;
    } else {
        q.mode = 1; q.s = s; q.r = 1.f / s;
    }
    return q;
}

// c = clamp(rne(w / s), qmin, qmax), decided on the exact quotient:
// k0 = rint(w * (1/s)) is within one of the answer; the signs of the exact
// residuals w - (k0 -+ 1/2) s (one fma each, exactly rounded, so the sign
// and zero-ness are exact) settle it, with ties to the even neighbour.
__device__ __forceinline__ int quant_code(float w, const QScale& q, int qmin, int qmax, int& bad) {
    if (q.mode == 0) { ++bad; return 0; }
    if (!(fabsf(w) <= 3.402823466e38f)) {
        ++bad;
        if (w != w) return 0;
        return w > 0.f ? qmax : qmin;
    }
    if (q.mode == 2) {
        if (fabsf(w) >= 0x1p60f) return w > 0.f ? qmax : qmin;  // |w/s| > 2^120
        w *= 0x1p64f;
    }
    float k0 = rintf(w * q.r);
    k0 = fminf(fmaxf(k0, (float)(qmin - 1)), (float)(qmax + 1));
    const float lo = fmaf(-(k0 - 0.5f), q.s, w);  // w - (k0 - 1/2) s
    const float hi = fmaf(-(k0 + 0.5f), q.s, w);  // w - (k0 + 1/2) s
    int k = (int)k0;
    const bool even = (k & 1) == 0;
    if (lo < 0.f) k -= 1;
    else if (lo == 0.f) k = even ? k : k - 1;
    else if (hi > 0.f) k += 1;
    else if (hi == 0.f) k = even ? k : k + 1;
    return min(max(k, qmin), qmax);
}

__device__ __forceinline__ void warp_count(int bad, int32_t* bad_count) {
    unsigned m = __activemask();
    int tot = bad;
#pragma unroll
    for (int o = 16; o; o >>= 1) tot += __shfl_xor_sync(m, tot, o);
    if (bad_count && (threadIdx.x & 31) == __ffs(m) - 1 && tot) atomicAdd(bad_count, tot);
}

// 2-bit container: one thread per uint32 word (16 codes).
template <int WT>
__global__ void __launch_bounds__(256) k_pack2(const void* __restrict__ W, int64_t N, int64_t K, int grid,
                                               const uint16_t* __restrict__ S, uint32_t* __restrict__ P,
                                               int32_t* __restrict__ bad_count) {
    const int64_t words_per_row = K / 16;
    const int64_t wi = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    int bad = 0;
    if (wi < N * words_per_row) {
        const int64_t n = wi / words_per_row, i = wi - n * words_per_row;
        const QScale q = make_qscale(S[n * (K / kGroup) + i / 8]);
        const int qmin = grid_qmin(grid), qmax = grid_qmax(grid), off = grid_offset(grid);
        uint32_t word = 0;
#pragma unroll
        for (int c4 = 0; c4 < 4; ++c4) {
            float v[4];
            WLoad<WT>::four(W, n * K + 16 * i + 4 * c4, v);
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const int k = 4 * c4 + e;  // code index in the word
                const uint32_t u = (uint32_t)(quant_code(v[e], q, qmin, qmax, bad) + off);
                word |= u << ((k & 1) ? 16 + (k - 1) : k);  // even -> bits 2m, odd -> bits 16+2m
            }
        }
        P[wi] = word;
    }
    warp_count(bad, bad_count);
}

// 3 bits: one thread per block of 32 codes (three bit-plane words).
template <int WT>
__global__ void __launch_bounds__(256) k_pack3(const void* __restrict__ W, int64_t N, int64_t K,
                                               const uint16_t* __restrict__ S, uint32_t* __restrict__ P,
                                               int32_t* __restrict__ bad_count) {
    const int64_t blocks_per_row = K / 32;
    const int64_t bi = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    int bad = 0;
    if (bi < N * blocks_per_row) {
        const int64_t n = bi / blocks_per_row, j = bi - n * blocks_per_row;
        const QScale q = make_qscale(S[n * (K / kGroup) + j / 4]);
        uint32_t p0 = 0, p1 = 0, p2 = 0;
#pragma unroll
        for (int c4 = 0; c4 < 8; ++c4) {
            float v[4];
            WLoad<WT>::four(W, n * K + 32 * j + 4 * c4, v);
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const int k = 4 * c4 + e;
                const uint32_t u = (uint32_t)(quant_code(v[e], q, -4, 3, bad) + 4);
                const int pos = (k & 1) ? 16 + (k >> 1) : (k >> 1);
                p0 |= (u & 1u) << pos;
                p1 |= ((u >> 1) & 1u) << pos;
                p2 |= ((u >> 2) & 1u) << pos;
            }
        }
        P[3 * bi + 0] = p0;
        P[3 * bi + 1] = p1;
        P[3 * bi + 2] = p2;
    }
    warp_count(bad, bad_count);
}

// 5 trits per byte (ternary): one thread per byte of the padded row.  Group
// byte b < 25 holds codes 5b .. 5b+4 of its group, byte 25 codes 125..127,
// as sum_i (c_i + 1) 3^i; padding bytes are written as zero.
template <int WT>
__global__ void __launch_bounds__(256) k_pack_b3(const void* __restrict__ W, int64_t N, int64_t K,
                                                 const uint16_t* __restrict__ S, uint8_t* __restrict__ P,
                                                 int32_t* __restrict__ bad_count) {
    const int64_t G = K / kGroup, RB = b3_row_bytes(K);
    const int64_t t = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    int bad = 0;
    if (t < N * RB) {
        const int64_t n = t / RB, a = t - n * RB;
        uint32_t v = 0;
        if (a < kB3GroupBytes * G) {
            const int64_t j = a / kB3GroupBytes;
            const int b = (int)(a - j * kB3GroupBytes);
            const QScale q = make_qscale(S[n * G + j]);
            const int64_t k0 = n * K + j * kGroup + 5 * b;
            uint32_t p3 = 1;
#pragma unroll
            for (int i = 0; i < 5; ++i) {
                if (i < 3 || b < 25) {
                    v += (uint32_t)(quant_code(WLoad<WT>::one(W, k0 + i), q, -1, 1, bad) + 1) * p3;
                    p3 *= 3u;
                }
            }
        }
        P[t] = (uint8_t)v;
    }
    warp_count(bad, bad_count);
}

// ---- unpack -------------------------------------------------------------------
__global__ void __launch_bounds__(256) k_unpack2(const uint32_t* __restrict__ P, int64_t nwords,
                                                 int8_t* __restrict__ C) {
    const int64_t wi = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (wi >= nwords) return;
    const uint32_t w = __ldg(P + wi);
    uint32_t out[4];
#pragma unroll
    for (int q = 0; q < 4; ++q) {
        uint32_t o = 0;
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            const int k = 4 * q + e;
            const int shift = (k & 1) ? 16 + (k - 1) : k;
            const int c = (int)((w >> shift) & 3u) - 2;
            o |= (uint32_t)(uint8_t)(int8_t)c << (8 * e);
        }
        out[q] = o;
    }
    reinterpret_cast<uint4*>(C)[wi] = make_uint4(out[0], out[1], out[2], out[3]);
}

__global__ void __launch_bounds__(256) k_unpack3(const uint32_t* __restrict__ P, int64_t nblocks,
                                                 int8_t* __restrict__ C) {
    const int64_t bi = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (bi >= nblocks) return;
    const uint32_t p0 = __ldg(P + 3 * bi), p1 = __ldg(P + 3 * bi + 1), p2 = __ldg(P + 3 * bi + 2);
    uint32_t out[8];
#pragma unroll
    for (int q = 0; q < 8; ++q) {
        uint32_t o = 0;
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            const int k = 4 * q + e;
            const int pos = (k & 1) ? 16 + (k >> 1) : (k >> 1);
            const uint32_t u = ((p0 >> pos) & 1u) | (((p1 >> pos) & 1u) << 1) | (((p2 >> pos) & 1u) << 2);
            o |= (uint32_t)(uint8_t)(int8_t)((int)u - 4) << (8 * e);
        }
        out[q] = o;
    }
    uint4* dst = reinterpret_cast<uint4*>(C) + 2 * bi;
    dst[0] = make_uint4(out[0], out[1], out[2], out[3]);
    dst[1] = make_uint4(out[4], out[5], out[6], out[7]);
}

// 5 trits per byte: one thread per group byte; digit i of byte value v is
// floor(v / 3^i) mod 3, the code that digit minus 1.
__global__ void __launch_bounds__(256) k_unpack_b3(const uint8_t* __restrict__ P, int64_t N, int64_t K,
                                                   int8_t* __restrict__ C) {
    const int64_t G = K / kGroup, RB = b3_row_bytes(K), per_row = kB3GroupBytes * G;
    const int64_t t = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (t >= N * per_row) return;
    const int64_t n = t / per_row, a = t - n * per_row;
    const int64_t j = a / kB3GroupBytes;
    const int b = (int)(a - j * kB3GroupBytes);
    uint32_t v = __ldg(P + n * RB + a);
    int8_t* out = C + n * K + j * kGroup + 5 * b;
#pragma unroll
    for (int i = 0; i < 5; ++i) {
        if (i < 3 || b < 25) {
            out[i] = (int8_t)((int)(v % 3u) - 1);
            v /= 3u;
        }
    }
}

inline unsigned nblk(int64_t threads) { return (unsigned)((threads + 255) / 256); }

}  // namespace

cudaError_t launch_scales(const void* W, int wt, int64_t N, int64_t K, int grid, uint16_t* S, cudaStream_t st) {
    const int64_t warps = N * (K / kGroup);
    const unsigned blocks = (unsigned)((warps + 7) / 8);
    if (wt == kF32) k_scales<kF32><<<blocks, 256, 0, st>>>(W, N, K, grid, S);
    else k_scales<kBF16><<<blocks, 256, 0, st>>>(W, N, K, grid, S);
    return cudaGetLastError();
}

cudaError_t launch_pack(const void* W, int wt, int64_t N, int64_t K, int grid, const uint16_t* S, void* P,
                        int32_t* bad_count, cudaStream_t st) {
    if (bad_count) {
        cudaError_t e = cudaMemsetAsync(bad_count, 0, sizeof(int32_t), st);
        if (e != cudaSuccess) return e;
    }
    uint32_t* out = static_cast<uint32_t*>(P);
    if (grid == kTernaryB3) {
        const int64_t n = N * b3_row_bytes(K);
        uint8_t* bytes = static_cast<uint8_t*>(P);
        if (wt == kF32) k_pack_b3<kF32><<<nblk(n), 256, 0, st>>>(W, N, K, S, bytes, bad_count);
        else k_pack_b3<kBF16><<<nblk(n), 256, 0, st>>>(W, N, K, S, bytes, bad_count);
    } else if (grid == kInt3) {
        const int64_t n = N * (K / 32);
        if (wt == kF32) k_pack3<kF32><<<nblk(n), 256, 0, st>>>(W, N, K, S, out, bad_count);
        else k_pack3<kBF16><<<nblk(n), 256, 0, st>>>(W, N, K, S, out, bad_count);
    } else {
        const int64_t n = N * (K / 16);
        if (wt == kF32) k_pack2<kF32><<<nblk(n), 256, 0, st>>>(W, N, K, grid, S, out, bad_count);
        else k_pack2<kBF16><<<nblk(n), 256, 0, st>>>(W, N, K, grid, S, out, bad_count);
    }
    return cudaGetLastError();
}

cudaError_t launch_unpack(const void* P, int grid, int64_t N, int64_t K, int8_t* C, cudaStream_t st) {
    const uint32_t* in = static_cast<const uint32_t*>(P);
    if (grid == kTernaryB3) {
        const int64_t n = N * kB3GroupBytes * (K / kGroup);
        k_unpack_b3<<<nblk(n), 256, 0, st>>>(static_cast<const uint8_t*>(P), N, K, C);
    } else if (grid == kInt3) {
        const int64_t n = N * (K / 32);
        k_unpack3<<<nblk(n), 256, 0, st>>>(in, n, C);
    } else {
        const int64_t n = N * (K / 16);
        k_unpack2<<<nblk(n), 256, 0, st>>>(in, n, C);
    }
    return cudaGetLastError();
}

}  // namespace tb
