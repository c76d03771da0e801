// tb_rowwarp.cu -- batch-1 GEMV in a single launch, one warp per output row:
// the 5-trits-per-byte ternary layout (every size), and the 2-bit container
// and 3-bit planes for problems small enough that the stream-K path's fixed
// cost (activation records, pipeline ramp, split-tile combine) would
// dominate.  y[n] = sum_j s[n][j] * sum_{k in group j} c[n][k] x[k].
//
// ThinkBit page "ThinkBit은 2비트 양자화에서 추론 능력 보존을 추론 평가로
// 검증한다" (onedev.kr/papers/1416), section 어떻게 동작하나: w = c * s, the
// per-layer grid, one bf16 scale per 128 weights.  The bit layouts are the
// library's (include/tb.h).
//
// One lane per 128-group (Z lanes per row, Z the smallest power of two >=
// the group count, at most 32; a warp serves 32 / Z rows at once when a row
// has fewer than 32 groups).  A lane reads its group's bytes (the warp's
// loads of one row are contiguous), turns each stored code u into the
// float c = u - offset exactly (2^23 + u as a float bit pattern, minus
// 2^23 + offset) and accumulates c * x in fp32 against the activations,
// which every CTA stages in shared memory as fp32, one padded row per
// group.  The group sum is scaled once; lanes of a row are combined by a
// fixed butterfly, so results are deterministic.
#include <algorithm>

#include "tb_device.cuh"
#include "tb_internal.h"

namespace tb {
namespace {

constexpr int kRWThreads = 256;
constexpr int kRWWarps = kRWThreads / 32;

// largest dynamic shared memory a CTA may use on sm_100a
constexpr size_t kRWMaxSmem = 227 * 1024;

// c = u - offset as a float, exact for small u
template <int OFF>
__device__ __forceinline__ float code_f(uint32_t u) {
    return __uint_as_float(0x4B000000u | u) - (8388608.0f + (float)OFF);
}

// One 128-group of one row: sum_k c_k x_k in fp32, k in order within each
// pair of codes the layout stores together.
template <int LAYOUT>
struct RowGroup;

// 5 trits per byte: 26 bytes, digit d = c + 1, byte b < 25 = codes 5b..5b+4,
// byte 25 = codes 125..127.  Staged rows of 129 floats: lanes on
// consecutive groups read consecutive banks with scalar loads.
template <>
struct RowGroup<kTernaryB3> {
    static constexpr int kStride = 129;
    static constexpr int kGroupBytes = (int)kB3GroupBytes;
    static __host__ __device__ int64_t row_bytes(int64_t K) { return b3_row_bytes(K); }
    static __device__ __forceinline__ float dot(const uint8_t* g, const float* xg) {
        // 26 j is even and rows start on 16 bytes: half-word loads are aligned
        const uint16_t* gp = reinterpret_cast<const uint16_t*>(g);
        float part = 0.f;
#pragma unroll
        for (int h = 0; h < 13; ++h) {
            const uint32_t w = __ldg(gp + h);  // group bytes 2h (low) and 2h + 1 (high)
#pragma unroll
            for (int e = 0; e < 2; ++e) {
                const int b = 2 * h + e;
                uint32_t v = e ? (w >> 8) : (w & 0xFFu);
#pragma unroll
                for (int i = 0; i < 5; ++i) {
                    if (i < 3 || b < 25) {                            // byte 25 holds three codes
                        const uint32_t q = __umulhi(v, 0x55555556u);  // floor(v / 3), v < 2^31
                        part = fmaf(code_f<1>(v - 3u * q), xg[5 * b + i], part);
                        v = q;
                    }
                }
            }
        }
        return part;
    }
};

// 2-bit container (ternary and 2-bit grids): 32 bytes = 8 words; in word q,
// code 16q+2m at bits 2m and code 16q+2m+1 at bits 16+2m: one shift and
// mask give both codes of the pair (k, k+1), read against x as a float2.
// Staged rows of 130 floats (8-byte aligned pairs; two wavefronts per load,
// the minimum for 64-bit loads).
template <>
struct RowGroup<kInt2> {
    static constexpr int kStride = 130;
    static constexpr int kGroupBytes = 32;
    static __host__ __device__ int64_t row_bytes(int64_t K) { return K / 4; }
    static __device__ __forceinline__ float dot(const uint8_t* g, const float* xg) {
        const uint4* p = reinterpret_cast<const uint4*>(g);  // 32 j: 16-byte aligned
        const uint4 a = __ldg(p), b = __ldg(p + 1);
        const uint32_t w[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
        float part = 0.f;
#pragma unroll
        for (int q = 0; q < 8; ++q) {
#pragma unroll
            for (int m = 0; m < 8; ++m) {
                const uint32_t t = (w[q] >> (2 * m)) & 0x00030003u;
                const float2 xv = *reinterpret_cast<const float2*>(xg + 16 * q + 2 * m);
                part = fmaf(code_f<2>(t & 0xFFFFu), xv.x, part);
                part = fmaf(code_f<2>(t >> 16), xv.y, part);
            }
        }
        return part;
    }
};

// 3 bits: 48 bytes = 4 blocks of planes p0 p1 p2; in block bq, code
// 32bq+2m is bit m of each plane and code 32bq+2m+1 bit 16+m.
template <>
struct RowGroup<kInt3> {
    static constexpr int kStride = 130;
    static constexpr int kGroupBytes = 48;
    static __host__ __device__ int64_t row_bytes(int64_t K) { return 3 * K / 8; }
    static __device__ __forceinline__ float dot(const uint8_t* g, const float* xg) {
        const uint4* p = reinterpret_cast<const uint4*>(g);  // 48 j: 16-byte aligned
        const uint4 a = __ldg(p), b = __ldg(p + 1), c = __ldg(p + 2);
        const uint32_t w[12] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w, c.x, c.y, c.z, c.w};
        float part = 0.f;
#pragma unroll
        for (int bq = 0; bq < 4; ++bq) {
            const uint32_t p0 = w[3 * bq], p1 = w[3 * bq + 1], p2 = w[3 * bq + 2];
#pragma unroll
            for (int m = 0; m < 16; ++m) {
                const uint32_t t = ((p0 >> m) & 0x00010001u) | (((p1 >> m) & 0x00010001u) << 1) |
                                   (((p2 >> m) & 0x00010001u) << 2);
                const float2 xv = *reinterpret_cast<const float2*>(xg + 32 * bq + 2 * m);
                part = fmaf(code_f<4>(t & 0xFFFFu), xv.x, part);
                part = fmaf(code_f<4>(t >> 16), xv.y, part);
            }
        }
        return part;
    }
};

template <int LAYOUT>
size_t rw_smem_bytes(int64_t K) {
    return (size_t)(K / kGroup) * RowGroup<LAYOUT>::kStride * sizeof(float);
}

template <int LAYOUT>
__global__ void __launch_bounds__(kRWThreads) k_gemv_rowwarp(const uint8_t* __restrict__ P,
                                                             const uint16_t* __restrict__ S,
                                                             const uint16_t* __restrict__ x, void* __restrict__ Y,
                                                             int ydt, int64_t N, int64_t K, int zlog) {
    constexpr int kStride = RowGroup<LAYOUT>::kStride;
    extern __shared__ __align__(16) float xs[];  // [G][kStride]
    const int G = (int)(K / kGroup);
    const int64_t RB = RowGroup<LAYOUT>::row_bytes(K);
    for (int64_t i = threadIdx.x; i < K; i += kRWThreads)
        xs[(i >> 7) * kStride + (i & 127)] = bf16_bits_to_float(__ldg(x + i));
    __syncthreads();

    const int lane = threadIdx.x & 31, Z = 1 << zlog, R = 32 >> zlog;
    const int r = lane >> zlog, jl = lane & (Z - 1);
    const int64_t wg = (int64_t)blockIdx.x * kRWWarps + (threadIdx.x >> 5);
    const int64_t stride = (int64_t)gridDim.x * kRWWarps * R;
    for (int64_t n0 = wg * R; n0 < N; n0 += stride) {  // warp-uniform
        const int64_t n = n0 + r;
        float acc = 0.f;
        if (n < N) {
            const uint8_t* row = P + n * RB;
            const uint16_t* srow = S + n * G;
            for (int j = jl; j < G; j += Z) {
                const float part = RowGroup<LAYOUT>::dot(row + RowGroup<LAYOUT>::kGroupBytes * j, xs + j * kStride);
                acc = fmaf(bf16_bits_to_float(__ldg(srow + j)), part, acc);
            }
        }
        for (int o = Z >> 1; o; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
        if (jl == 0 && n < N) {
            if (ydt == kF32) static_cast<float*>(Y)[n] = acc;
            else static_cast<__nv_bfloat16*>(Y)[n] = __float2bfloat16_rn(acc);
        }
    }
}

template <int LAYOUT>
cudaError_t launch_rowwarp(const void* packed, const uint16_t* scales, const uint16_t* x, void* y, int ydt, int64_t N,
                           int64_t K, cudaStream_t st) {
    static bool ready[64] = {false};
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
    if (!ready[dev]) {
        e = cudaFuncSetAttribute((const void*)k_gemv_rowwarp<LAYOUT>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 (int)kRWMaxSmem);
        if (e != cudaSuccess) return e;
        ready[dev] = true;
    }
    const size_t smem = rw_smem_bytes<LAYOUT>(K);
    const int64_t G = K / kGroup;
    int zlog = 0;
    while ((1 << zlog) < G && zlog < 5) ++zlog;
    const int64_t rows_per_warp_step = 32 >> zlog;
    int sms = 0, per_sm = 0;
    if ((e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess) return e;
    if ((e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, k_gemv_rowwarp<LAYOUT>, kRWThreads, smem)) !=
        cudaSuccess)
        return e;
    if (per_sm < 1) return cudaErrorInvalidConfiguration;
    const int64_t want = (N + kRWWarps * rows_per_warp_step - 1) / (kRWWarps * rows_per_warp_step);
    const int64_t ctas = std::max<int64_t>(1, std::min<int64_t>(want, (int64_t)sms * per_sm));
    k_gemv_rowwarp<LAYOUT><<<(unsigned)ctas, kRWThreads, smem, st>>>(static_cast<const uint8_t*>(packed), scales, x,
                                                                       y, ydt, N, K, zlog);
    return cudaGetLastError();
}

}  // namespace

bool gemv_rowwarp_supported(int grid, int64_t K) {
    switch (grid) {
        case kTernaryB3: return rw_smem_bytes<kTernaryB3>(K) <= kRWMaxSmem;
        case kInt3: return rw_smem_bytes<kInt3>(K) <= kRWMaxSmem;
        default: return rw_smem_bytes<kInt2>(K) <= kRWMaxSmem;
    }
}

cudaError_t launch_gemv_rowwarp(const void* packed, int grid, const uint16_t* scales, const uint16_t* x, void* y,
                                int ydt, int64_t N, int64_t K, cudaStream_t st) {
    switch (grid) {
        case kTernaryB3: return launch_rowwarp<kTernaryB3>(packed, scales, x, y, ydt, N, K, st);
        case kInt3: return launch_rowwarp<kInt3>(packed, scales, x, y, ydt, N, K, st);
        default: return launch_rowwarp<kInt2>(packed, scales, x, y, ydt, N, K, st);  // ternary and 2-bit
    }
}

}  // namespace tb
